"""Pins of the CPU oracle against what the pages and the mathematics fix.

Each pin is chosen so that a plausible slip in the oracle (a dropped term, a
wrong sign, group or centroid index, a transposed operand, a wrong bit order)
fails at least one test:

* packing: hand-derived golden rows (bit order, nibble order, 3-bit word
  straddles) and round trips;
* Eq. 1 (SpaLLM, section 2.2): fancy-index dequantisation equals the literal
  one-hot sketching matrix product, and Pi has exactly one 1 per row;
* the identity example (SpaLLM, section 2.4): a full-rank identity held
  exactly by the two shared values {0, 1};
* a dense special case (group size = k, idx[i, j] = j mod k) that reduces every
  product to a library matmul;
* the corrected Eq. 6 ("Sketch to Adapt" discussion, reply Q1): the binned
  gradient equals dY (M X)^T computed through M, obeys the partition
  invariant, and equals central finite differences of L = sum(Y * dY);
* task routing (SpaLLM, section 2.3): LUT sets are independent per token;
* the counts the pages print (22M trainables, 160M LoRA, >= 32x).
"""
import os

import numpy as np
import pytest

import oracle
from compressive_fine_tuning_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# ---------------------------------------------------------------------------
# packing
# ---------------------------------------------------------------------------

def _read_pack_fixtures():
    rows = []
    with open(os.path.join(GOLDEN, "pack_layout.txt")) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            bits, d, spec, hexbytes = [p.strip() for p in line.split("|")]
            bits, d = int(bits), int(d)
            idx = np.zeros(d, dtype=np.uint8)
            if spec == "ramp16":
                idx[:] = np.arange(d) % 16
            elif spec == "ramp4":
                idx[:] = np.arange(d) % 4
            else:
                for item in spec.split():
                    j, v = item.split(":")
                    idx[int(j)] = int(v)
            expect = np.array([int(h, 16) for h in hexbytes.split()], dtype=np.uint8)
            rows.append((bits, d, idx, expect))
    return rows


PACK_FIXTURES = _read_pack_fixtures()


@pytest.mark.parametrize("bits,d,idx,expect", PACK_FIXTURES)
def test_pack_golden(bits, d, idx, expect):
    got = oracle.pack(idx[None, :], bits)
    assert got.shape == (1, expect.size)
    np.testing.assert_array_equal(got[0], expect)
    np.testing.assert_array_equal(oracle.unpack(expect[None, :], 1, d, bits)[0], idx)


def test_pack_fixture_count():
    assert len(PACK_FIXTURES) == 5
    assert {b for b, *_ in PACK_FIXTURES} == {2, 3, 4}


@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("d", [32, 96, 160, 1376])
def test_pack_roundtrip(bits, d):
    rng = synth.rng_for(100 + bits + d)
    idx = rng.integers(0, 1 << bits, size=(5, d), dtype=np.uint8)
    p = oracle.pack(idx, bits)
    assert p.shape == (5, oracle.row_stride_bytes(d, bits))
    assert p.shape[1] % 16 == 0
    np.testing.assert_array_equal(oracle.unpack(p, 5, d, bits), idx)
    # the padding past the data is zero
    used = (d * bits + 7) // 8
    assert not p[:, used:].any()


def test_pack_every_3bit_straddle():
    # each index alone at its maximum value, one row per position
    idx = np.zeros((32, 64), dtype=np.uint8)
    for j in range(32):
        idx[j, j] = 7
        idx[j, 32 + (31 - j)] = 5
    p = oracle.pack(idx, 3)
    np.testing.assert_array_equal(oracle.unpack(p, 32, 64, 3), idx)
    # three set bits per lone 7, two per lone 5
    assert all(int(np.unpackbits(p[j]).sum()) == 5 for j in range(32))


def test_row_stride():
    assert oracle.row_stride_bytes(4096, 4) == 2048
    assert oracle.row_stride_bytes(11008, 4) == 5504
    assert oracle.row_stride_bytes(11008, 2) == 2752
    assert oracle.row_stride_bytes(5120, 3) == 1920
    assert oracle.row_stride_bytes(13824, 3) == 5184
    assert oracle.row_stride_bytes(96, 2) == 32      # 24 data bytes padded to 32
    assert oracle.row_stride_bytes(32, 3) == 16      # 12 data bytes padded to 16


# ---------------------------------------------------------------------------
# Eq. 1 with groups per row
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("gpr", [1, 2, 4])
@pytest.mark.parametrize("bits", [2, 3, 4])
def test_dequant_is_pi_times_w(gpr, bits):
    c = synth.layer_case(7, n=6, d=64, bits=bits, gpr=gpr, T=1)
    a = oracle.dequant(c.idx, c.lut[0])
    b = oracle.dequant_via_sketch_matrix(c.idx, c.lut[0])
    np.testing.assert_array_equal(a, b)


def test_sketch_matrix_one_hot_rows():
    c = synth.layer_case(8, n=4, d=64, bits=4, gpr=2, T=1)
    gs = 32
    for i in range(4):
        for g in range(2):
            pi = oracle.sketch_matrix(c.idx[i, g * gs:(g + 1) * gs], 16)
            assert pi.shape == (gs, 16)
            np.testing.assert_array_equal(pi.sum(axis=1), np.ones(gs))
            assert set(np.unique(pi)) <= {0.0, 1.0}
    cnt = oracle.bin_counts(c.idx, 2, 16)
    np.testing.assert_array_equal(cnt.sum(axis=2), np.full((4, 2), gs))


def test_dequant_group_boundary():
    # columns 0..15 use group 0's table and 16..31 group 1's, nothing else
    idx = np.zeros((1, 32), dtype=np.uint8)
    lut = np.zeros((1, 2, 4), dtype=np.float16)
    lut[0, 0, 0] = 1.0
    lut[0, 1, 0] = -2.0
    th = oracle.dequant(idx, lut)
    np.testing.assert_array_equal(th[0, :16], 1.0)
    np.testing.assert_array_equal(th[0, 16:], -2.0)


# ---------------------------------------------------------------------------
# identity example (SpaLLM, section 2.4)
# ---------------------------------------------------------------------------

def identity_case(n, T, seed=3):
    rng = synth.rng_for(seed)
    idx = np.eye(n, dtype=np.uint8)            # 1 on the diagonal, 0 elsewhere
    lut = np.full((1, n, 1, 4), np.nan, dtype=np.float16)
    lut[..., 0] = 0.0
    lut[..., 1] = 1.0                            # entries 2, 3 are never selected
    x = synth.bf16_bits_to_f64(synth.make_bf16(rng, (T, n), 1.0))
    dy = synth.bf16_bits_to_f64(synth.make_bf16(rng, (T, n), 1e-2))
    return idx, lut, x, dy


@pytest.mark.parametrize("n", [64, 512])
def test_identity_two_values(n):
    idx, lut, x, dy = identity_case(n, T=5)
    np.testing.assert_array_equal(oracle.dequant(idx, lut[0]), np.eye(n))
    np.testing.assert_array_equal(oracle.forward(x, idx, lut), x)
    np.testing.assert_array_equal(oracle.backward_input(dy, idx, lut), dy)
    dw = oracle.backward_lut(x, dy, idx, 1, 4)
    np.testing.assert_allclose(dw[:, 0, 1], (dy * x).sum(axis=0), rtol=1e-12, atol=0)
    total = dy.T @ x
    np.testing.assert_allclose(dw[:, 0, 0], total.sum(axis=1) - np.diag(total), rtol=1e-9, atol=1e-12)
    np.testing.assert_array_equal(dw[:, 0, 2:], 0.0)


# ---------------------------------------------------------------------------
# dense special case: group size = k and idx[i, j] = j mod k lays the LUT out
# as an arbitrary dense matrix, so every product is a library matmul
# ---------------------------------------------------------------------------

def dense_case(n=24, d=64, T=7, ntask=1, seed=11):
    rng = synth.rng_for(seed)
    k = 16
    gpr = d // k
    idx = np.tile(np.arange(d) % k, (n, 1)).astype(np.uint8)
    lut = rng.normal(0, 0.05, size=(ntask, n, gpr, k)).astype(np.float16)
    x = synth.bf16_bits_to_f64(synth.make_bf16(rng, (T, d), 1.0))
    dy = synth.bf16_bits_to_f64(synth.make_bf16(rng, (T, n), 1e-2))
    return idx, lut, x, dy, gpr, k


def test_dense_forward_is_matmul():
    idx, lut, x, dy, gpr, k = dense_case()
    theta = lut[0].astype(np.float64).reshape(idx.shape)   # [n, d]
    np.testing.assert_allclose(oracle.forward(x, idx, lut), np.matmul(x, theta.T), rtol=1e-12, atol=1e-14)


def test_dense_backward_input_is_matmul():
    idx, lut, x, dy, gpr, k = dense_case()
    theta = lut[0].astype(np.float64).reshape(idx.shape)
    np.testing.assert_allclose(oracle.backward_input(dy, idx, lut), np.matmul(dy, theta), rtol=1e-12, atol=1e-16)


def test_dense_backward_lut_is_dense_gradient():
    idx, lut, x, dy, gpr, k = dense_case()
    dw = oracle.backward_lut(x, dy, idx, gpr, k)
    np.testing.assert_allclose(dw.reshape(idx.shape), np.matmul(dy.T, x), rtol=1e-12, atol=1e-16)


# ---------------------------------------------------------------------------
# the corrected Eq. 6
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("gpr,bits", [(1, 2), (2, 3), (4, 4)])
def test_eq6_routes_agree(gpr, bits):
    c = synth.layer_case(21, n=10, d=64, bits=bits, gpr=gpr, T=6)
    np.testing.assert_allclose(oracle.eq6_forward(c.x, c.idx, c.lut[0]),
                               oracle.forward(c.x, c.idx, c.lut), rtol=1e-12, atol=1e-15)
    np.testing.assert_allclose(oracle.eq6_backward_lut(c.x, c.dy, c.idx, gpr, c.k),
                               oracle.backward_lut(c.x, c.dy, c.idx, gpr, c.k), rtol=1e-10, atol=1e-15)


@pytest.mark.parametrize("gpr", [1, 2])
def test_partition_invariant(gpr):
    c = synth.layer_case(22, n=12, d=128, bits=3, gpr=gpr, T=9)
    dw = oracle.backward_lut(c.x, c.dy, c.idx, gpr, c.k)
    dense = np.matmul(c.dy.T, c.x).reshape(12, gpr, 128 // gpr).sum(axis=2)
    np.testing.assert_allclose(dw.sum(axis=2), dense, rtol=1e-10, atol=1e-14)


def _loss(x, idx, lut, dy, task=None):
    return float((oracle.forward(x, idx, lut, task) * dy).sum())


def test_lut_gradient_finite_differences():
    c = synth.layer_case(23, n=5, d=64, bits=2, gpr=2, T=4)
    lut = c.lut.astype(np.float64)
    dw = oracle.backward_lut(c.x, c.dy, c.idx, c.gpr, c.k)
    h = 1e-3
    fd = np.zeros_like(dw)
    for i in range(c.n):
        for g in range(c.gpr):
            for cc in range(c.k):
                lp = lut.copy(); lp[0, i, g, cc] += h
                lm = lut.copy(); lm[0, i, g, cc] -= h
                fd[i, g, cc] = (_loss(c.x, c.idx, lp, c.dy) - _loss(c.x, c.idx, lm, c.dy)) / (2 * h)
    # L is linear in w, so central differences are exact up to rounding
    np.testing.assert_allclose(fd, dw, rtol=1e-7, atol=1e-11)


def test_input_gradient_finite_differences():
    c = synth.layer_case(24, n=6, d=32, bits=4, gpr=1, T=3)
    dx = oracle.backward_input(c.dy, c.idx, c.lut)
    h = 1e-3
    fd = np.zeros_like(dx)
    for t in range(c.T):
        for j in range(c.d):
            xp = c.x.copy(); xp[t, j] += h
            xm = c.x.copy(); xm[t, j] -= h
            fd[t, j] = (_loss(xp, c.idx, c.lut, c.dy) - _loss(xm, c.idx, c.lut, c.dy)) / (2 * h)
    np.testing.assert_allclose(fd, dx, rtol=1e-7, atol=1e-12)


def test_lut_gradient_sign_and_scale():
    # one token, one row, one column: dw[0, 0, idx] = dy * x exactly
    idx = np.array([[2] + [0] * 31], dtype=np.uint8)
    x = np.zeros((1, 32)); x[0, 0] = 3.0
    dy = np.array([[-0.5]])
    dw = oracle.backward_lut(x, dy, idx, 1, 4)
    expect = np.zeros((1, 1, 4)); expect[0, 0, 2] = -1.5
    np.testing.assert_array_equal(dw, expect)


# ---------------------------------------------------------------------------
# several LUT sets sharing one index map (SpaLLM, section 2.3)
# ---------------------------------------------------------------------------

def test_task_routing_is_per_token():
    c = synth.layer_case(31, n=8, d=64, bits=4, gpr=2, T=10, ntask=3)
    y = oracle.forward(c.x, c.idx, c.lut, c.task)
    dx = oracle.backward_input(c.dy, c.idx, c.lut, c.task)
    for t in range(c.T):
        tau = int(c.task[t])
        one = c.lut[tau:tau + 1]
        np.testing.assert_allclose(y[t], oracle.forward(c.x[t:t + 1], c.idx, one)[0], rtol=1e-13, atol=0)
        np.testing.assert_allclose(dx[t], oracle.backward_input(c.dy[t:t + 1], c.idx, one)[0], rtol=1e-13, atol=0)
    dw = oracle.backward_lut(c.x, c.dy, c.idx, c.gpr, c.k, task=c.task, ntask=3)
    for tau in range(3):
        rows = c.task == tau
        np.testing.assert_allclose(dw[tau], oracle.backward_lut(c.x[rows], c.dy[rows], c.idx, c.gpr, c.k),
                                   rtol=1e-12, atol=1e-15)


def test_task_ids_validated():
    c = synth.layer_case(32, n=4, d=32, bits=2, gpr=1, T=3, ntask=2)
    with pytest.raises(ValueError):
        oracle.forward(c.x, c.idx, c.lut, np.array([0, 2, 1], dtype=np.int32))
    with pytest.raises(ValueError):
        oracle.forward(c.x, c.idx, c.lut, None)


# ---------------------------------------------------------------------------
# counts printed on the pages
# ---------------------------------------------------------------------------

def _read_counts():
    out = {}
    with open(os.path.join(GOLDEN, "paper_counts.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                p = [s.strip() for s in line.split("|")]
                out[p[0]] = (float(p[5]), float(p[6]))
    return out


def test_page_counts():
    counts = _read_counts()
    v, tol = counts["spallm_gpr1_4bit_trainables"]
    got = oracle.trainable_params(synth.LLAMA2_7B, 32, 1, 16)
    assert got == 21_757_952 and abs(got - v) <= tol
    v, tol = counts["lora_r64_trainables"]
    got = oracle.lora_params(synth.LLAMA2_7B, 32, 64)
    assert got == 159_907_840 and abs(got - v) <= tol
    v, _ = counts["min_compression_factor_7b"]
    factors = [oracle.compression_factor(c, g, k) for c in (4096, 11008) for g in (1, 2, 4, 8) for k in (4, 8, 16)]
    assert min(factors) == v
    v, tol = counts["llama3_70b_4bit_gpr4_bytes"]
    got = oracle.sketched_model_bytes(synth.LLAMA3_70B, 80, 4, 4, dense_params=2 * 128256 * 8192)
    idx_bytes = 80 * sum(n * d for n, d in synth.LLAMA3_70B) // 2
    assert idx_bytes == 34_225_520_640 and abs(got - v) <= tol


# ---------------------------------------------------------------------------
# the input recipe itself
# ---------------------------------------------------------------------------

def test_synth_recipe():
    for bits in (2, 3, 4):
        b = synth.base_lut(bits).astype(np.float64)
        assert b.size == 1 << bits and np.all(np.diff(b) > 0)
        np.testing.assert_allclose(b, -b[::-1], rtol=0, atol=0)   # symmetric quantiles
    cent = np.array([-1.0, 0.0, 2.0], dtype=np.float16)
    got = synth.nearest_centroid(np.array([-0.5, -0.4, 1.0, 1.01, 5.0, -9.0]), cent)
    np.testing.assert_array_equal(got, [0, 1, 1, 2, 2, 0])          # ties go low
    bits16 = synth.f32_to_bf16_bits(np.array([1.0, 1.00390625, 1.01171875, -2.0], dtype=np.float32))
    np.testing.assert_array_equal(bits16, [0x3F80, 0x3F80, 0x3F82, 0xC000])  # RNE
