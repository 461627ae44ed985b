"""Helpers shared by the GPU parity tests: move seeded cases to the device,
and the tolerance checks (fp32 accumulation, bf16 weights and bf16 outputs)."""
from __future__ import annotations

import numpy as np
import torch

import oracle
from compressive_fine_tuning_b200 import synth

# Y and dX: the per-element bound  |err| <= 1e-2 * ||ref row||_2  and a tighter
# gate  |err| <= 2^-8 * (|X| |Theta_hat|^T) + 2^-8 * |ref|  that covers the bf16
# rounding of each weight (relative 2^-9) and of the output (2^-9) with a
# factor-two margin; fp32 accumulation error is orders of magnitude smaller.
ROW_TOL = 1e-2
GATE = 2.0 ** -8
# dlut: ||err||_F <= 2e-3 ||ref||_F and, per (row, group),
# ||err||_2 <= 2e-3 ||ref[i, g]||_2 + 1e-6 ||ref||_inf
DLUT_REL = 2e-3


def dev_case(c: synth.LayerCase, device="cuda"):
    from compressive_fine_tuning_b200 import sk
    idx = torch.from_numpy(c.idx).to(device)
    packed = sk.pack(idx, c.bits)
    lut = torch.from_numpy(c.lut).to(device)
    X = torch.from_numpy(c.x_bits.view(np.int16)).to(device).view(torch.bfloat16)
    dY = torch.from_numpy(c.dy_bits.view(np.int16)).to(device).view(torch.bfloat16)
    task = None if c.task is None else torch.from_numpy(c.task).to(device)
    return packed, lut, X, dY, task


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    bits = t.detach().contiguous().view(torch.int16).cpu().numpy().view(np.uint16)
    return synth.bf16_bits_to_f64(bits)


def check_rows(got: np.ndarray, ref: np.ndarray, absbound: np.ndarray, what: str):
    err = np.abs(got - ref)
    row = np.linalg.norm(ref, axis=1, keepdims=True)
    bad = err > ROW_TOL * row + 1e-30
    assert not bad.any(), f"{what}: {bad.sum()} elements beyond 1e-2*||row||; worst {err.max():.3e}"
    gate = GATE * absbound + GATE * np.abs(ref) + 1e-30
    bad = err > gate
    assert not bad.any(), (f"{what}: {bad.sum()} elements beyond the bf16 gate; "
                           f"worst ratio {(err / gate).max():.3f} at {np.unravel_index((err / gate).argmax(), err.shape)}")


def check_fwd(c: synth.LayerCase, Y: torch.Tensor, rows=None):
    idx, lut = c.idx, c.lut
    if rows is not None:
        idx, lut = idx[rows], lut[:, rows]
    ref = oracle.forward(c.x, idx, lut, c.task)
    bound = oracle.forward(np.abs(c.x), idx, np.abs(lut.astype(np.float64)), c.task)
    got = bf16_to_f64(Y)
    if rows is not None:
        got = got[:, rows]
    check_rows(got, ref, bound, "Y")


def check_bwd_input(c: synth.LayerCase, dX: torch.Tensor):
    ref = oracle.backward_input(c.dy, c.idx, c.lut, c.task)
    bound = oracle.backward_input(np.abs(c.dy), c.idx, np.abs(c.lut.astype(np.float64)), c.task)
    check_rows(bf16_to_f64(dX), ref, bound, "dX")


def check_dlut(got: np.ndarray, ref: np.ndarray, what="dlut"):
    got = np.asarray(got, dtype=np.float64).reshape(ref.shape)
    fro = np.linalg.norm(ref)
    err = np.linalg.norm(got - ref)
    assert err <= DLUT_REL * fro + 1e-30, f"{what}: relative Frobenius error {err / max(fro, 1e-300):.3e}"
    per = np.linalg.norm(got - ref, axis=-1)
    lim = DLUT_REL * np.linalg.norm(ref, axis=-1) + 1e-6 * np.abs(ref).max()
    bad = per > lim
    assert not bad.any(), f"{what}: {bad.sum()} (row, group) bins beyond tolerance"
