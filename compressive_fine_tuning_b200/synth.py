"""Seeded synthetic inputs for the sketched linear layer.

This module only draws inputs.  It holds none of the layer's arithmetic (no
dequantisation, no matmul, no binning), so both the CPU oracle under
``oracle/`` and the CUDA path can be fed from it without sharing any of the
method.

Recipe (restating the workloads of "SpaLLM: Unified Compressive Adaptation of
LLMs with Sketching", section 2.2 and section 3, on LLaMA-shaped layers):

* base LUT: the ``k = 2**bits`` centroids are sorted Gaussian quantiles
  ``0.02 * Phi^-1((c + 0.5) / k)``, computed in float64 and rounded to fp16
  (round-to-nearest-even);
* index map: ``theta ~ N(0, 0.02)`` drawn in float64 and mapped to the nearest
  base centroid (ties to the lowest centroid), which stands in for the
  sketching stage that the pages run on real weights;
* per-(task, row, group) LUTs: the base LUT times a seeded factor
  ``U(0.5, 1.5)`` rounded to fp16, a stand-in for fine-tuned tables (identical
  tables would hide row, group and task indexing mistakes);
* activations ``X ~ N(0, 1)`` and output gradients ``dY ~ N(0, 0.01)``
  (second parameter = standard deviation), rounded to bf16;
* task ids uniform over ``[0, ntask)``.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np
from scipy.special import ndtri

LUT_STD = 0.02
X_STD = 1.0
DY_STD = 1e-2


def rng_for(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round-to-nearest-even); return raw uint16 bits."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    u = x.view(np.uint32)
    # u + 0x7FFF + (bit 16 of u), in uint32: finite inputs stay below 2^32
    # (the largest finite pattern is 0xFF7FFFFF)
    t = u >> np.uint32(16)
    t &= np.uint32(1)
    t += np.uint32(0x7FFF)
    t += u
    t >>= np.uint32(16)
    r = t.astype(np.uint16)
    nan = np.isnan(x)
    if nan.any():
        r[nan] = 0x7FC0
    return r


def bf16_bits_to_f64(b: np.ndarray) -> np.ndarray:
    """Widen raw bf16 bits exactly to float64."""
    u = (np.asarray(b, dtype=np.uint16).astype(np.uint32) << 16)
    return u.view(np.float32).astype(np.float64)


def base_lut(bits: int, std: float = LUT_STD) -> np.ndarray:
    """Sorted Gaussian-quantile centroids, fp16, shape [k]."""
    k = 1 << bits
    q = ndtri((np.arange(k, dtype=np.float64) + 0.5) / k) * std
    return q.astype(np.float16)


def nearest_centroid(theta: np.ndarray, centroids_f16: np.ndarray) -> np.ndarray:
    """Index of the nearest centroid for each theta (ties to the lowest index).

    ``centroids_f16`` must be sorted ascending and distinct.  A value exactly on
    a midpoint goes to the lower centroid: the answer is the number of
    midpoints strictly below theta.
    """
    v = centroids_f16.astype(np.float64)
    assert np.all(np.diff(v) > 0)
    mid = (v[:-1] + v[1:]) * 0.5  # exact in float64 for fp16 inputs
    return np.searchsorted(mid, theta, side="left").astype(np.uint8)


def make_idx(rng: np.random.Generator, n: int, d: int, bits: int,
             chunk_rows: int = 1024) -> np.ndarray:
    """uint8 [n, d] index map: nearest base centroid of theta ~ N(0, 0.02)."""
    cent = base_lut(bits)
    out = np.empty((n, d), dtype=np.uint8)
    for r0 in range(0, n, chunk_rows):
        r1 = min(n, r0 + chunk_rows)
        theta = rng.normal(0.0, LUT_STD, size=(r1 - r0, d))
        out[r0:r1] = nearest_centroid(theta, cent)
    return out


def make_lut(rng: np.random.Generator, ntask: int, n: int, gpr: int, bits: int,
             jitter: bool = True) -> np.ndarray:
    """fp16 [ntask, n, gpr, k] LUTs: base centroids times a seeded U(0.5, 1.5) factor."""
    base = base_lut(bits).astype(np.float64)
    if not jitter:
        return np.broadcast_to(base.astype(np.float16), (ntask, n, gpr, base.size)).copy()
    f = rng.uniform(0.5, 1.5, size=(ntask, n, gpr, 1))
    return (f * base[None, None, None, :]).astype(np.float16)


def make_bf16(rng: np.random.Generator, shape, std: float) -> np.ndarray:
    """Raw bf16 bits (uint16) of N(0, std) samples."""
    return f32_to_bf16_bits(rng.normal(0.0, std, size=shape).astype(np.float32))


def make_task(rng: np.random.Generator, T: int, ntask: int) -> np.ndarray:
    return rng.integers(0, ntask, size=T, dtype=np.int32)


@dataclasses.dataclass
class LayerCase:
    """One sketched linear layer and one batch of activations / gradients."""
    n: int
    d: int
    bits: int
    gpr: int
    T: int
    ntask: int
    idx: np.ndarray            # uint8 [n, d]
    lut: np.ndarray            # fp16 [ntask, n, gpr, k]
    x_bits: np.ndarray         # uint16 (bf16) [T, d]
    dy_bits: np.ndarray        # uint16 (bf16) [T, n]
    task: Optional[np.ndarray]  # int32 [T] or None (single LUT set)

    @property
    def k(self) -> int:
        return 1 << self.bits

    @property
    def x(self) -> np.ndarray:
        return bf16_bits_to_f64(self.x_bits)

    @property
    def dy(self) -> np.ndarray:
        return bf16_bits_to_f64(self.dy_bits)


def layer_case(seed: int, n: int, d: int, bits: int, gpr: int, T: int,
               ntask: int = 1, jitter: bool = True, with_task: Optional[bool] = None) -> LayerCase:
    rng = rng_for(seed)
    idx = make_idx(rng, n, d, bits)
    lut = make_lut(rng, ntask, n, gpr, bits, jitter=jitter)
    x = make_bf16(rng, (T, d), X_STD)
    dy = make_bf16(rng, (T, n), DY_STD)
    if with_task is None:
        with_task = ntask > 1
    task = make_task(rng, T, ntask) if with_task else None
    return LayerCase(n, d, bits, gpr, T, ntask, idx, lut, x, dy, task)


# LLaMA-shaped layer lists (n = out features, d = in features).
LLAMA2_7B = [(4096, 4096)] * 4 + [(11008, 4096)] * 2 + [(4096, 11008)]
LLAMA2_13B = [(5120, 5120)] * 4 + [(13824, 5120)] * 2 + [(5120, 13824)]
LLAMA3_70B = [(8192, 8192), (1024, 8192), (1024, 8192), (8192, 8192),
              (28672, 8192), (28672, 8192), (8192, 28672)]
LAYER_NAMES = ["q_proj", "k_proj", "v_proj", "o_proj", "gate_proj", "up_proj", "down_proj"]


# ---------------------------------------------------------------------------
# Sketching-stage inputs ("SpaLLM", section 2.2: dense weights and a small
# calibration set of layer inputs; the pages use 128 sequences of 2048 tokens)
# ---------------------------------------------------------------------------

CALIB_COL_SIGMA = 0.5


@dataclasses.dataclass
class SketchCase:
    """A dense weight and calibration activations for the sketching stage."""
    n: int
    d: int
    s: int
    theta: np.ndarray       # float32 [n, d], N(0, 0.02)
    x_bits: np.ndarray      # uint16 (bf16) [s, d]

    @property
    def x(self) -> np.ndarray:
        return bf16_bits_to_f64(self.x_bits)


def make_calib(rng: np.random.Generator, s: int, d: int) -> np.ndarray:
    """Raw bf16 bits [s, d]: N(0, 1) activations times a per-column scale
    exp(N(0, 0.5)), so that columns differ in energy as layer inputs do."""
    scale = np.exp(rng.normal(0.0, CALIB_COL_SIGMA, size=(1, d)))
    return f32_to_bf16_bits((rng.normal(0.0, 1.0, size=(s, d)) * scale).astype(np.float32))


def sketch_case(seed: int, n: int, d: int, s: int) -> SketchCase:
    rng = rng_for(seed)
    theta = rng.normal(0.0, LUT_STD, size=(n, d)).astype(np.float32)
    return SketchCase(n, d, s, theta, make_calib(rng, s, d))


def make_upper(rng: np.random.Generator, d: int) -> np.ndarray:
    """float64 [d, d] upper-triangular matrix with a positive diagonal
    (U(0.5, 1.5)) and N(0, 0.3 / sqrt(d)) entries above it: an arbitrary
    inverse-Hessian factor for testing the mapping step on its own."""
    u = np.triu(rng.normal(0.0, 0.3 / np.sqrt(d), size=(d, d)), 1)
    u[np.diag_indices(d)] = rng.uniform(0.5, 1.5, size=d)
    return u


def make_hinv_diag(rng: np.random.Generator, d: int) -> np.ndarray:
    """float64 [d] positive inverse-Hessian diagonals spread over two decades."""
    return 10.0 ** rng.uniform(-1.0, 1.0, size=d)
