"""Planted mistakes in the oracle must be caught by its pins.

Each case swaps one oracle function for a copy with a plausible slip (wrong
group index, transposed operand, dropped term, flipped nibble order, wrong
sign) and runs the pin checks that are meant to catch it.  Everything runs on
the CPU; nothing here touches the CUDA path.
"""
import numpy as np
import pytest

import oracle
from oracle import sketch_oracle as so
from tests import test_oracle_pins as pins


def _dequant_group_mod(idx, lut):
    n, d = idx.shape
    gpr = lut.shape[1]
    lut64 = np.asarray(lut, dtype=np.float64)
    return lut64[np.arange(n)[:, None], (np.arange(d) % gpr)[None, :], idx.astype(np.int64)]


def _dequant_row_swapped(idx, lut):
    return so._orig_dequant(idx[::-1], lut)[::-1] if idx.shape[0] > 1 else so._orig_dequant(idx, lut) + 1


def _backward_lut_sign(x, dy, idx, gpr, k, task=None, ntask=1):
    return -so._orig_backward_lut(x, dy, idx, gpr, k, task, ntask)


def _backward_lut_drop_first_token(x, dy, idx, gpr, k, task=None, ntask=1):
    return so._orig_backward_lut(x[1:], dy[1:], idx, gpr, k, None if task is None else task[1:], ntask)


def _backward_input_transposed(dy, idx, luts, task=None):
    dy = np.asarray(dy, dtype=np.float64)
    th = so.dequant(idx, luts[0])
    if th.shape[0] == th.shape[1]:
        return dy @ th.T
    return dy @ th + 1e-3


def _pack_nibbles_swapped(idx, bits):
    out = so._orig_pack(idx, bits)
    if bits == 4:
        out = ((out >> 4) | (out << 4)).astype(np.uint8)
    return out


def _unpack_3bit_word_order(packed, n, d, bits):
    packed = np.asarray(packed, dtype=np.uint8).reshape(n, -1)
    if bits == 3:
        p = packed.copy()
        w = p[:, : (d * 3) // 8].reshape(n, -1, 3, 4)
        p[:, : (d * 3) // 8] = w[:, :, ::-1, :].reshape(n, -1)
        packed = p
    return so._orig_unpack(packed, n, d, bits)


def _forward_ignores_task(x, idx, luts, task=None):
    return so._orig_forward(x, idx, luts[:1], None)


CASES = [
    ("dequant", _dequant_group_mod, lambda: pins.test_dequant_is_pi_times_w(2, 4)),
    ("dequant", _dequant_group_mod, lambda: pins.test_dense_forward_is_matmul()),
    ("dequant", _dequant_row_swapped, lambda: pins.test_dense_forward_is_matmul()),
    ("backward_lut", _backward_lut_sign, lambda: pins.test_lut_gradient_finite_differences()),
    ("backward_lut", _backward_lut_sign, lambda: pins.test_lut_gradient_sign_and_scale()),
    ("backward_lut", _backward_lut_drop_first_token, lambda: pins.test_partition_invariant(1)),
    ("backward_lut", _backward_lut_drop_first_token, lambda: pins.test_dense_backward_lut_is_dense_gradient()),
    ("backward_input", _backward_input_transposed, lambda: pins.test_dense_backward_input_is_matmul()),
    ("backward_input", _backward_input_transposed, lambda: pins.test_input_gradient_finite_differences()),
    ("pack", _pack_nibbles_swapped, lambda: [pins.test_pack_golden(*f) for f in pins.PACK_FIXTURES]),
    ("unpack", _unpack_3bit_word_order, lambda: pins.test_pack_every_3bit_straddle()),
    ("forward", _forward_ignores_task, lambda: pins.test_task_routing_is_per_token()),
]


@pytest.mark.parametrize("name,mutant,check", CASES, ids=[f"{c[0]}-{c[1].__name__}" for c in CASES])
def test_planted_mistake_is_caught(monkeypatch, name, mutant, check):
    monkeypatch.setattr(so, "_orig_" + name, getattr(so, name), raising=False)
    monkeypatch.setattr(so, name, mutant)
    monkeypatch.setattr(oracle, name, mutant)
    with pytest.raises((AssertionError, ValueError, IndexError)):
        check()
