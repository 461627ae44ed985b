"""Parity of the LUT update kernels (bin counts, AdamW, SGD) with the oracle.

Bin counts are integers and must match bit for bit.  The updates run in fp32
on the device and in fp64 in the oracle: master values and moments must agree
to a few fp32 ulps over several steps, and the fp16 LUTs the layer reads to
within one fp16 ulp (the fp32 master may sit on the other side of an fp16
rounding tie).
"""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

import oracle  # noqa: E402
from compressive_fine_tuning_b200 import synth  # noqa: E402
from tests import gpu_cases as gc  # noqa: E402

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from compressive_fine_tuning_b200 import sk  # noqa: F401
    yield
    torch.cuda.synchronize()


@pytest.mark.parametrize("bits,n,d,gpr", [(2, 8, 64, 1), (3, 40, 1376, 43), (4, 136, 320, 5), (4, 64, 4096, 8)])
def test_bin_counts_exact(bits, n, d, gpr):
    from compressive_fine_tuning_b200 import sk
    c = synth.layer_case(42000 + bits + n, n=n, d=d, bits=bits, gpr=gpr, T=1)
    packed, *_ = gc.dev_case(c)
    got = sk.bin_counts(packed, bits, gpr, n, d).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.bin_counts(c.idx, gpr, 1 << bits))
    assert (got.sum(axis=-1) == d // gpr).all()


def _close(got, want, what):
    np.testing.assert_allclose(got, want, rtol=2e-5, atol=1e-6 * (np.abs(want).max() + 1e-30), err_msg=what)


def _fp16_within_one_ulp(lut16, master64):
    """Every fp16 LUT value is within one fp16 spacing of the oracle's value."""
    a = np.asarray(lut16, dtype=np.float16).astype(np.float64)
    b = np.asarray(master64, dtype=np.float64).astype(np.float16).astype(np.float64)
    tol = np.spacing(np.maximum(np.abs(a), np.abs(b)).astype(np.float16)).astype(np.float64)
    assert (np.abs(a - b) <= tol).all(), float(np.max(np.abs(a - b) - tol))


@pytest.mark.parametrize("averaged", [False, True])
@pytest.mark.parametrize("wd", [0.0, 0.01])
def test_adamw_matches_oracle(averaged, wd):
    from compressive_fine_tuning_b200 import sk
    bits, ntask, n, d, gpr = 4, 2, 48, 512, 4
    c = synth.layer_case(42100, n=n, d=d, bits=bits, gpr=gpr, T=1)
    packed, *_ = gc.dev_case(c)
    counts = sk.bin_counts(packed, bits, gpr, n, d) if averaged else None
    counts_np = oracle.bin_counts(c.idx, gpr, 16) if averaged else None
    rng = synth.rng_for(42101)
    shape = (ntask, n, gpr, 16)
    p = (rng.standard_normal(shape) * 0.02 + 0.2).astype(np.float32)
    master = torch.from_numpy(p.copy()).cuda()
    m = torch.zeros_like(master)
    v = torch.zeros_like(master)
    lut = torch.empty(shape, dtype=torch.float16, device="cuda")
    P, M, V = p.astype(np.float64), np.zeros(shape), np.zeros(shape)
    lr, b1, b2, eps = 1e-3, 0.9, 0.99, 1e-8
    for step in range(1, 4):
        g = (rng.standard_normal(shape) * 1e-3).astype(np.float32)
        sk.lut_adamw_(master, m, v, torch.from_numpy(g).cuda(), bits, step, lr, b1, b2, eps, wd, counts=counts, lut=lut)
        P, M, V = oracle.adamw_step(P, M, V, g, step, lr, b1, b2, eps, wd, counts=counts_np)
        _close(master.cpu().numpy(), P, "master")
        _close(m.cpu().numpy(), M, "m")
        _close(v.cpu().numpy(), V, "v")
        _fp16_within_one_ulp(lut.cpu().numpy(), P)


def test_sgd_matches_oracle():
    from compressive_fine_tuning_b200 import sk
    bits, n, gpr = 2, 16, 2
    rng = synth.rng_for(42200)
    shape = (3, n, gpr, 4)
    p = (rng.standard_normal(shape) * 0.1).astype(np.float32)
    g = (rng.standard_normal(shape)).astype(np.float32)
    master = torch.from_numpy(p.copy()).cuda()
    lut = torch.empty(shape, dtype=torch.float16, device="cuda")
    sk.lut_sgd_(master, torch.from_numpy(g).cuda(), bits, 0.01, lut=lut)
    want = oracle.sgd_step(p, g, 0.01)
    _close(master.cpu().numpy(), want, "master")
    _fp16_within_one_ulp(lut.cpu().numpy(), want)


def test_one_training_step_end_to_end():
    """forward -> loss sum(Y * dY) -> LUT gradient -> AdamW -> forward again,
    on the device and in the oracle; the second forward must meet the usual
    Y bounds against the oracle's updated LUTs."""
    from compressive_fine_tuning_b200 import sk
    c = synth.layer_case(42300, n=256, d=1024, bits=4, gpr=4, T=96)
    packed, lut16, X, dY, task = gc.dev_case(c)
    master = lut16.float().contiguous()
    m, v = torch.zeros_like(master), torch.zeros_like(master)
    grad = sk.linear_bwd_lut(packed, 4, 4, X, dY, None, 1)
    sk.lut_adamw_(master, m, v, grad.reshape(master.shape).contiguous(), 4, 1, 1e-3, lut=lut16)
    # oracle: the same step in fp64 from the same fp16 LUT, then rounded to fp16
    g_ref = oracle.backward_lut(c.x, c.dy, c.idx, 4, 16)[None]
    P, _, _ = oracle.adamw_step(c.lut.astype(np.float64), np.zeros(g_ref.shape), np.zeros(g_ref.shape), g_ref, 1,
                                1e-3, 0.9, 0.999, 1e-8, 0.0)
    new_lut = lut16.cpu().numpy()
    _fp16_within_one_ulp(new_lut, P)
    c2 = synth.LayerCase(c.n, c.d, c.bits, c.gpr, c.T, c.ntask, c.idx, new_lut, c.x_bits, c.dy_bits, None)
    gc.check_fwd(c2, sk.linear_fwd(packed, lut16, 4, X, None))
