"""Parity of the sketching-stage kernels with the oracle (SpaLLM section 2.2).

* Gram matrix: fp32 tensor-core accumulation of s products against the
  float64 oracle, per element within s * 2^-23 * sqrt(H_ii H_jj): the
  worst-case bound of fp32 summation (unit roundoff 2^-23 covers an
  accumulator that truncates) times sum_t |x_ti x_tj| <= sqrt(H_ii H_jj).
* Inverse factor: float64 on both sides from the same fp32 H; U and
  diag(H^-1) within 1e-9 relative to their largest entries.
* Lloyd and the mapping make integer decisions against float32 midpoints and
  carry float64 sums on both sides, so LUTs (fp16 bits), update counts and
  index maps must match exactly given the same inputs.
* The whole chain with the GPU's own Gram matrix differs from the oracle's
  float64 Gram matrix in the last fp32 bits, so it is checked by properties:
  almost all LUT entries and indices identical, and the same output error.
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from compressive_fine_tuning_b200 import synth  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from compressive_fine_tuning_b200 import sk  # noqa: F401
    yield
    torch.cuda.synchronize()


def _sk():
    from compressive_fine_tuning_b200 import sk
    return sk


def _bf16(bits_u16: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(bits_u16.view(np.int16)).cuda().view(torch.bfloat16)


def _check_word():
    return _sk().device_check(clear=True)


# ---------------------------------------------------------------------------
# Gram matrix
# ---------------------------------------------------------------------------

def _check_gram(got: np.ndarray, want: np.ndarray, s: int):
    dg = np.sqrt(np.abs(np.diag(want)))
    bound = s * 2.0 ** -23 * dg[:, None] * dg[None, :] + 1e-30
    err = np.abs(got - want)
    assert (err <= bound).all(), f"worst ratio {(err / bound).max():.3f}"


@pytest.mark.parametrize("s,d", [(1, 64), (64, 64), (1000, 136), (777, 520), (4100, 1024)])
def test_gram_matches_oracle(s, d):
    c = synth.make_calib(synth.rng_for(60000 + s + d), s, d)
    H = _sk().gram(_bf16(c))
    _check_gram(H.cpu().double().numpy(), oracle.gram(synth.bf16_bits_to_f64(c)), s)
    assert _check_word() == 0


def test_gram_accumulates_batches():
    rng = synth.rng_for(60001)
    a, b = synth.make_calib(rng, 300, 192), synth.make_calib(rng, 517, 192)
    H = _sk().gram(_bf16(a))
    _sk().gram(_bf16(b), H, accumulate=True)
    want = oracle.gram(synth.bf16_bits_to_f64(np.concatenate([a, b])))
    _check_gram(H.cpu().double().numpy(), want, 817)


def test_gram_of_no_tokens():
    X = torch.empty((0, 128), dtype=torch.bfloat16, device="cuda")
    H = torch.full((128, 128), 7.0, device="cuda")
    _sk().gram(X, H, accumulate=True)
    assert (H == 7.0).all()
    _sk().gram(X, H)
    assert (H == 0.0).all()


def test_gram_full_size_sampled():
    """The calibration set of the pages (128 x 2048 tokens) on a 4096-wide
    layer input; 96 sampled entries against float64 dot products."""
    s, d = 128 * 2048, 4096
    g = torch.Generator(device="cuda").manual_seed(60002)
    X = torch.randn((s, d), generator=g, device="cuda", dtype=torch.float32).to(torch.bfloat16)
    H = _sk().gram(X)
    rng = synth.rng_for(60003)
    ii, jj = rng.integers(0, d, 96), rng.integers(0, d, 96)
    ii[:8] = jj[:8]                                           # a few diagonal entries
    Xi = X[:, torch.from_numpy(ii).cuda()].double()
    Xj = X[:, torch.from_numpy(jj).cuda()].double()
    want = (Xi * Xj).sum(0).cpu().numpy()
    got = H[torch.from_numpy(ii).cuda(), torch.from_numpy(jj).cuda()].double().cpu().numpy()
    dg = X.float().pow(2).sum(0).double().cpu().numpy()
    bound = s * 2.0 ** -23 * np.sqrt(dg[ii] * dg[jj])
    assert (np.abs(got - want) <= bound).all()
    del X, H
    torch.cuda.empty_cache()


# ---------------------------------------------------------------------------
# Inverse factor
# ---------------------------------------------------------------------------

def _gram_f32(seed, d, s=None):
    x = synth.bf16_bits_to_f64(synth.make_calib(synth.rng_for(seed), s or 3 * d, d))
    return oracle.gram(x).astype(np.float32)


@pytest.mark.parametrize("d", [1, 40, 64, 65, 200, 331, 1024])
def test_inverse_factor_matches_oracle(d):
    h32 = _gram_f32(60010 + d, d)
    U, hd = _sk().inverse_factor(torch.from_numpy(h32).cuda(), 0.01)
    u_ref, hd_ref = oracle.inverse_factor(oracle.damped(np.triu(h32.astype(np.float64)) +
                                                        np.triu(h32.astype(np.float64), 1).T, 0.01))
    U = U.cpu().numpy()
    assert np.all(np.tril(U, -1) == 0.0)
    np.testing.assert_allclose(U, u_ref, rtol=0, atol=1e-9 * np.abs(u_ref).max())
    np.testing.assert_allclose(hd.cpu().numpy(), hd_ref, rtol=1e-9)
    assert _check_word() == 0


def test_inverse_factor_dead_column_and_upper_triangle_only():
    d = 96
    h = _gram_f32(60020, d).astype(np.float64)
    h[:, 17] = 0.0
    h[17, :] = 0.0
    h_in = np.triu(h) + np.tril(np.full((d, d), np.nan), -1)    # the lower triangle is never read
    U, hd = _sk().inverse_factor(torch.from_numpy(h_in.astype(np.float32)).cuda(), 0.05)
    u_ref, hd_ref = oracle.inverse_factor(oracle.damped(h, 0.05))
    np.testing.assert_allclose(U.cpu().numpy(), u_ref, rtol=0, atol=1e-9 * np.abs(u_ref).max())
    np.testing.assert_allclose(hd.cpu().numpy(), hd_ref, rtol=1e-9)


def test_inverse_factor_flags_a_matrix_that_is_not_positive_definite():
    h = -np.eye(64, dtype=np.float32)
    _sk().inverse_factor(torch.from_numpy(h).cuda(), 0.0)
    assert _check_word() & _sk().SK_CHECK_NOT_SPD


def test_inverse_factor_full_size():
    """A 4096-wide layer input: the factor of the damped fp32 Gram matrix."""
    d = 4096
    h32 = _gram_f32(60030, d, 2 * d)
    U, hd = _sk().inverse_factor(torch.from_numpy(h32).cuda(), 0.01)
    h = h32.astype(np.float64)
    u_ref, hd_ref = oracle.inverse_factor(oracle.damped(np.triu(h) + np.triu(h, 1).T, 0.01))
    np.testing.assert_allclose(U.cpu().numpy(), u_ref, rtol=0, atol=1e-8 * np.abs(u_ref).max())
    np.testing.assert_allclose(hd.cpu().numpy(), hd_ref, rtol=1e-8)
    assert _check_word() == 0


# ---------------------------------------------------------------------------
# Weighted Lloyd
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits,n,d,gpr", [(2, 8, 64, 1), (3, 12, 96, 1), (4, 24, 1024, 8), (4, 10, 1376, 1),
                                          (2, 6, 4096, 2), (3, 3, 2000, 5)])
def test_lloyd_matches_oracle(bits, n, d, gpr):
    rng = synth.rng_for(60100 + bits * 7 + d)
    theta = (rng.standard_normal((n, d)) * 0.02).astype(np.float32)
    hd = synth.make_hinv_diag(rng, d)
    lut, iters = _sk().lloyd(torch.from_numpy(theta).cuda(), torch.from_numpy(hd).cuda(), bits, gpr, 100)
    want = oracle.lloyd_luts(theta, hd, bits, gpr, 100)
    np.testing.assert_array_equal(lut.cpu().numpy().view(np.uint16), want.view(np.uint16))
    gs = d // gpr
    it_ref = [[oracle.lloyd(theta[i, g * gs:(g + 1) * gs], hd[g * gs:(g + 1) * gs], 1 << bits, 100)[2]
               for g in range(gpr)] for i in range(n)]
    np.testing.assert_array_equal(iters.cpu().numpy(), np.array(it_ref))


@pytest.mark.parametrize("max_iter", [0, 1, 3])
def test_lloyd_iteration_cap(max_iter):
    rng = synth.rng_for(60200 + max_iter)
    theta = (rng.standard_normal((5, 512)) * 0.02).astype(np.float32)
    hd = synth.make_hinv_diag(rng, 512)
    lut, iters = _sk().lloyd(torch.from_numpy(theta).cuda(), torch.from_numpy(hd).cuda(), 4, 2, max_iter)
    want = oracle.lloyd_luts(theta, hd, 4, 2, max_iter)
    np.testing.assert_array_equal(lut.cpu().numpy().view(np.uint16), want.view(np.uint16))
    assert (iters.cpu().numpy() <= max_iter).all()


def test_lloyd_longest_group_and_constant_groups():
    rng = synth.rng_for(60300)
    theta = (rng.standard_normal((3, 16384)) * 0.02).astype(np.float32)
    theta[2] = 0.0125                                  # a constant row
    hd = synth.make_hinv_diag(rng, 16384)
    lut, _ = _sk().lloyd(torch.from_numpy(theta).cuda(), torch.from_numpy(hd).cuda(), 4, 1, 100)
    want = oracle.lloyd_luts(theta, hd, 4, 1, 100)
    np.testing.assert_array_equal(lut.cpu().numpy().view(np.uint16), want.view(np.uint16))


def test_lloyd_full_size_sampled():
    """Every group of a 4096 x 4096 layer (GPR = 8, 4-bit); 48 sampled groups
    against the oracle."""
    n, d, gpr, bits = 4096, 4096, 8, 4
    rng = synth.rng_for(60400)
    theta = (rng.standard_normal((n, d)) * 0.02).astype(np.float32)
    hd = synth.make_hinv_diag(rng, d)
    lut, iters = _sk().lloyd(torch.from_numpy(theta).cuda(), torch.from_numpy(hd).cuda(), bits, gpr, 100)
    lut = lut.cpu().numpy().view(np.uint16)
    gs = d // gpr
    for e in rng.integers(0, n * gpr, 48):
        i, g = divmod(int(e), gpr)
        cent, _, _ = oracle.lloyd(theta[i, g * gs:(g + 1) * gs], hd[g * gs:(g + 1) * gs], 1 << bits, 100)
        np.testing.assert_array_equal(lut[i, g], cent.astype(np.float16).view(np.uint16))


# ---------------------------------------------------------------------------
# Mapping with error compensation
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits,n,d,gpr", [(2, 5, 32, 1), (4, 40, 200, 5), (3, 17, 256, 2), (4, 64, 1024, 8),
                                          (2, 33, 520, 4), (3, 7, 195, 3), (4, 129, 65, 1)])
def test_sketch_round_matches_oracle(bits, n, d, gpr):
    rng = synth.rng_for(60500 + n + d)
    theta = (rng.standard_normal((n, d)) * 0.02).astype(np.float32)
    u = synth.make_upper(rng, d)
    lut = synth.make_lut(rng, 1, n, gpr, bits)[0]
    idx = _sk().sketch_round(torch.from_numpy(theta).cuda(), torch.from_numpy(u).cuda(),
                             torch.from_numpy(lut).cuda(), bits)
    np.testing.assert_array_equal(idx.cpu().numpy(), oracle.sketch_round(theta, u, lut))
    assert _check_word() == 0


def test_sketch_round_flags_a_descending_lut():
    rng = synth.rng_for(60600)
    theta = (rng.standard_normal((4, 64)) * 0.02).astype(np.float32)
    lut = synth.make_lut(rng, 1, 4, 1, 2)[0][..., ::-1].copy()
    _sk().sketch_round(torch.from_numpy(theta).cuda(), torch.from_numpy(np.eye(64)).cuda(),
                       torch.from_numpy(lut).cuda(), 2)
    assert _check_word() & _sk().SK_CHECK_LUT_ORDER


def test_sketch_round_full_size_sampled_rows():
    """A 4096 x 4096 layer; rows are independent given U and their LUTs, so
    16 sampled rows are mapped by the oracle and compared."""
    n, d, gpr, bits = 4096, 4096, 8, 4
    rng = synth.rng_for(60700)
    theta = (rng.standard_normal((n, d)) * 0.02).astype(np.float32)
    u = synth.make_upper(rng, d)
    lut = synth.make_lut(rng, 1, n, gpr, bits)[0]
    idx = _sk().sketch_round(torch.from_numpy(theta).cuda(), torch.from_numpy(u).cuda(),
                             torch.from_numpy(lut).cuda(), bits).cpu().numpy()
    rows = rng.choice(n, 16, replace=False)
    np.testing.assert_array_equal(idx[rows], oracle.sketch_round(theta[rows], u, lut[rows]))


# ---------------------------------------------------------------------------
# The whole stage
# ---------------------------------------------------------------------------

def test_chain_from_a_shared_gram_matrix_matches_exactly():
    """inverse factor -> Lloyd -> mapping on the device from the same fp32 H
    the oracle uses: LUTs and index map identical."""
    n, d, gpr, bits = 48, 512, 4, 4
    c = synth.sketch_case(60800, n, d, 2048)
    h32 = oracle.gram(c.x).astype(np.float32)
    packed, lut, idx = _sk().sketch_layer(torch.from_numpy(c.theta).cuda(), None, bits, gpr,
                                          H=torch.from_numpy(h32).cuda())
    u_ref, hd_ref = oracle.inverse_factor(oracle.damped(h32.astype(np.float64), 0.01))
    lut_ref = oracle.lloyd_luts(c.theta, hd_ref, bits, gpr, 100)
    idx_ref = oracle.sketch_round(c.theta, u_ref, lut_ref)
    np.testing.assert_array_equal(lut.cpu().numpy().view(np.uint16), lut_ref.view(np.uint16))
    np.testing.assert_array_equal(idx.cpu().numpy(), idx_ref)
    np.testing.assert_array_equal(packed.cpu().numpy(), oracle.pack(idx_ref, bits))


def test_chain_with_device_gram_matches_by_properties():
    n, d, gpr, bits = 64, 512, 2, 3
    c = synth.sketch_case(60900, n, d, 4096)
    _, lut, idx = _sk().sketch_layer(torch.from_numpy(c.theta).cuda(), _bf16(c.x_bits), bits, gpr)
    idx_ref, lut_ref = oracle.sketch_layer(c.theta, c.x, bits, gpr)
    lut, idx = lut.cpu().numpy(), idx.cpu().numpy()
    assert (lut == lut_ref).mean() >= 0.99
    assert (idx == idx_ref).mean() >= 0.98
    h = oracle.damped(oracle.gram(c.x), 0.01)
    got = oracle.proxy_loss(c.theta, oracle.dequant(idx, lut), h)
    want = oracle.proxy_loss(c.theta, oracle.dequant(idx_ref, lut_ref), h)
    assert abs(got - want) <= 0.01 * want


@pytest.mark.parametrize("bits", [2, 4])
def test_identity_is_sketched_exactly_on_the_device(bits):
    """SpaLLM section 2.4: the identity is represented exactly by two values."""
    d = 128
    x = synth.make_calib(synth.rng_for(61000), 512, d)
    packed, lut, idx = _sk().sketch_layer(torch.eye(d, device="cuda"), _bf16(x), bits, 1)
    np.testing.assert_array_equal(oracle.dequant(idx.cpu().numpy(), lut.cpu().numpy()), np.eye(d))


def test_sketched_linear_module_from_dense():
    """SketchedLinear.from_dense runs the stage on the device; its forward and
    LUT gradient match the oracle evaluated on the module's own index map and
    LUTs, two LUT sets route per token, and the gradient of the fp32 master
    LUTs is the unrounded fp32 LUT gradient (dY ~ N(0, 1e-2), 1024 tokens,
    the 2e-3 bounds of the parity tests)."""
    from tests import gpu_cases as gc
    sk = _sk()
    n, d, gpr, bits, T = 128, 256, 2, 4, 1024
    c = synth.sketch_case(61100, n, d, 1024)
    mod = sk.SketchedLinear.from_dense(torch.from_numpy(c.theta).cuda(), _bf16(c.x_bits), bits, gpr, ntask=2)
    assert mod.lut.dtype == torch.float32 and mod.lut16.dtype == torch.float16
    idx = sk.unpack(mod.packed, n, d, bits).cpu().numpy()
    lut = mod.lut16.cpu().numpy()
    np.testing.assert_array_equal(mod.lut.detach().cpu().numpy(), lut.astype(np.float32))
    rng = synth.rng_for(61101)
    xb = synth.make_bf16(rng, (T, d), synth.X_STD)
    dyb = synth.make_bf16(rng, (T, n), synth.DY_STD)
    task = synth.make_task(rng, T, 2)
    X = _bf16(xb)
    Y = mod(X, torch.from_numpy(task).cuda())
    x64 = synth.bf16_bits_to_f64(xb)
    ref = oracle.forward(x64, idx, lut, task)
    absb = oracle.forward(np.abs(x64), idx, np.abs(lut.astype(np.float64)), task)
    gc.check_rows(gc.bf16_to_f64(Y), ref, absb, "module forward")
    Y.backward(_bf16(dyb))
    assert mod.lut.grad.dtype == torch.float32
    dl_ref = oracle.backward_lut(x64, synth.bf16_bits_to_f64(dyb), idx, gpr, 1 << bits, task=task, ntask=2)
    gc.check_dlut(mod.lut.grad.cpu().numpy(), dl_ref, "module lut.grad (fp32)")

    # a torch optimizer changes the master in place: the fp16 tables follow it
    with torch.no_grad():
        mod.lut.mul_(1.25)
    Y2 = mod(X, torch.from_numpy(task).cuda())
    lut2 = mod.lut16.cpu().numpy()
    np.testing.assert_array_equal(lut2, (mod.lut.detach().cpu().numpy()).astype(np.float16))
    gc.check_rows(gc.bf16_to_f64(Y2), oracle.forward(x64, idx, lut2, task),
                  oracle.forward(np.abs(x64), idx, np.abs(lut2.astype(np.float64)), task), "module forward after step")
    # the library's AdamW step rewrites master and fp16 tables together
    m, v = torch.zeros_like(mod.lut), torch.zeros_like(mod.lut)
    mod.adamw_step(m, v, step=1, lr=1e-3)
    np.testing.assert_array_equal(mod.lut16.cpu().numpy(), mod.lut.detach().cpu().numpy().astype(np.float16))
