"""Parity of the CUDA path (through the C ABI) with the CPU oracle.

Integer work (pack, unpack, dequantised bf16 weights) must match bit for bit;
Y and dX must meet the per-row bound and the bf16 gate in gpu_cases; the LUT
gradient must meet the 2e-3 relative bounds.  Shapes span several tiles with
ragged tails; token counts cross every dispatch threshold.
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
    from compressive_fine_tuning_b200 import sk  # noqa: F401  (fails loudly if the library is missing)
    torch.manual_seed(0)
    yield
    torch.cuda.synchronize()


def _sk():
    from compressive_fine_tuning_b200 import sk
    return sk


# ---------------------------------------------------------------------------
# a0 / a1: packing and dequantisation, bit-exact
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 3, 4])
@pytest.mark.parametrize("n,d", [(1, 32), (37, 96), (40, 1376), (9, 4096)])
def test_pack_unpack_bit_exact(bits, n, d):
    sk = _sk()
    rng = synth.rng_for(1000 + 7 * bits + d)
    idx = rng.integers(0, 1 << bits, size=(n, d), dtype=np.uint8)
    got = sk.pack(torch.from_numpy(idx).cuda(), bits).cpu().numpy()
    np.testing.assert_array_equal(got, oracle.pack(idx, bits))
    back = sk.unpack(torch.from_numpy(oracle.pack(idx, bits)).cuda(), n, d, bits).cpu().numpy()
    np.testing.assert_array_equal(back, idx)
    assert sk.device_check() == 0


def test_pack_flags_out_of_range_index():
    sk = _sk()
    idx = np.zeros((8, 64), dtype=np.uint8)
    idx[3, 5] = 17   # 4-bit index out of range
    sk.device_check(clear=True)
    got = sk.pack(torch.from_numpy(idx).cuda(), 4).cpu().numpy()
    assert sk.device_check(clear=True) & sk.SK_CHECK_INDEX_RANGE
    masked = idx.copy(); masked[3, 5] = 17 & 15
    np.testing.assert_array_equal(got, oracle.pack(masked, 4))


@pytest.mark.parametrize("bits,gpr", [(2, 1), (2, 8), (3, 1), (3, 4), (4, 1), (4, 8), (4, 43)])
def test_dequant_bit_exact(bits, gpr):
    sk = _sk()
    d = 1376 if gpr == 43 else 512
    if gpr == 8 and d % (32 * gpr):
        d = 2048
    c = synth.layer_case(2000 + bits * 10 + gpr, n=48, d=d, bits=bits, gpr=gpr, T=1, ntask=2)
    packed, lut, *_ = gc.dev_case(c)
    for task in (0, 1):
        got = sk.dequant(packed, lut, bits, c.d, task).view(torch.int16).cpu().numpy().view(np.uint16)
        ref = synth.f32_to_bf16_bits(oracle.dequant(c.idx, c.lut[task]).astype(np.float32))
        np.testing.assert_array_equal(got, ref)


# ---------------------------------------------------------------------------
# a2-a4: forward, input gradient, LUT gradient
# ---------------------------------------------------------------------------

SHAPES = [
    # n, d, bits, gpr
    (256, 512, 4, 1),      # the tiny configuration
    (136, 320, 2, 5),      # ragged n and d, 64-column groups
    (264, 1376, 3, 1),     # one 1376-column group (down_proj-like group size)
    (128, 2752, 4, 2),     # 1376-column groups, two per row
    (64, 512, 4, 16),      # 32-column groups
    (200, 640, 2, 2),
]
TOKENS = [1, 3, 16, 67, 300]


def _case(shape, T, seed, ntask=1):
    n, d, bits, gpr = shape
    return synth.layer_case(seed, n=n, d=d, bits=bits, gpr=gpr, T=T, ntask=ntask)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("T", TOKENS)
def test_forward(shape, T):
    sk = _sk()
    c = _case(shape, T, 3000 + T)
    packed, lut, X, dY, task = gc.dev_case(c)
    Y = sk.linear_fwd(packed, lut, c.bits, X, task)
    gc.check_fwd(c, Y)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("T", TOKENS)
def test_bwd_input(shape, T):
    sk = _sk()
    c = _case(shape, T, 4000 + T)
    packed, lut, X, dY, task = gc.dev_case(c)
    dX = sk.linear_bwd_input(packed, lut, c.bits, c.d, dY, task)
    gc.check_bwd_input(c, dX)


@pytest.mark.parametrize("shape", SHAPES)
@pytest.mark.parametrize("T", TOKENS)
def test_bwd_lut(shape, T):
    sk = _sk()
    c = _case(shape, T, 5000 + T)
    packed, lut, X, dY, task = gc.dev_case(c)
    dl = sk.linear_bwd_lut(packed, c.bits, c.gpr, X, dY, task, 1)
    ref = oracle.backward_lut(c.x, c.dy, c.idx, c.gpr, c.k)
    gc.check_dlut(dl.cpu().numpy()[0], ref)


def test_bwd_lut_accumulate():
    sk = _sk()
    c = _case((128, 512, 4, 2), 20, 5100)
    packed, lut, X, dY, task = gc.dev_case(c)
    base = torch.full((1, c.n, c.gpr, c.k), 0.25, dtype=torch.float32, device="cuda")
    sk.linear_bwd_lut(packed, c.bits, c.gpr, X, dY, None, 1, out=base, accumulate=True)
    ref = oracle.backward_lut(c.x, c.dy, c.idx, c.gpr, c.k) + 0.25
    gc.check_dlut(base.cpu().numpy()[0], ref)


# ---------------------------------------------------------------------------
# several LUT sets (SpaLLM section 2.3)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("T", [1, 7, 64, 300])
def test_multitask(T):
    sk = _sk()
    c = synth.layer_case(6000 + T, n=128, d=1024, bits=4, gpr=4, T=T, ntask=8)
    packed, lut, X, dY, task = gc.dev_case(c)
    gc.check_fwd(c, sk.linear_fwd(packed, lut, c.bits, X, task))
    gc.check_bwd_input(c, sk.linear_bwd_input(packed, lut, c.bits, c.d, dY, task))
    dl = sk.linear_bwd_lut(packed, c.bits, c.gpr, X, dY, task, 8)
    ref = oracle.backward_lut(c.x, c.dy, c.idx, c.gpr, c.k, task=c.task, ntask=8)
    gc.check_dlut(dl.cpu().numpy(), ref)
    assert sk.device_check() == 0


def test_task_id_out_of_range_is_flagged():
    sk = _sk()
    c = synth.layer_case(6100, n=64, d=256, bits=4, gpr=1, T=5, ntask=3)
    c.task[2] = 7
    packed, lut, X, dY, task = gc.dev_case(c)
    sk.device_check(clear=True)
    Y = sk.linear_fwd(packed, lut, c.bits, X, task)
    assert sk.device_check(clear=True) & sk.SK_CHECK_TASK_RANGE
    assert float(Y[2].abs().max()) == 0.0
    ok = np.array([0, 1, 3, 4])
    sub = synth.LayerCase(c.n, c.d, c.bits, c.gpr, 4, c.ntask, c.idx, c.lut, c.x_bits[ok], c.dy_bits[ok], c.task[ok])
    gc.check_fwd(sub, Y[torch.from_numpy(ok).cuda()])


# ---------------------------------------------------------------------------
# pinned special cases
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n", [512, 4096])
@pytest.mark.parametrize("T", [1, 16, 300])
def test_identity_exact(n, T):
    """SpaLLM section 2.4: the identity held by two shared values is exact,
    so Y == X and dX == dY bit for bit (the unused entries are NaN)."""
    sk = _sk()
    rng = synth.rng_for(7000 + n + T)
    idx = torch.eye(n, dtype=torch.uint8, device="cuda")
    packed = sk.pack(idx, 2)
    lut = torch.full((1, n, 1, 4), float("nan"), dtype=torch.float16, device="cuda")
    lut[..., 0] = 0.0
    lut[..., 1] = 1.0
    X = torch.from_numpy(synth.make_bf16(rng, (T, n), 1.0).view(np.int16)).cuda().view(torch.bfloat16)
    dY = torch.from_numpy(synth.make_bf16(rng, (T, n), 1e-2).view(np.int16)).cuda().view(torch.bfloat16)
    Y = sk.linear_fwd(packed, lut, 2, X)
    assert torch.equal(Y.view(torch.int16), X.view(torch.int16))
    dX = sk.linear_bwd_input(packed, lut, 2, n, dY)
    assert torch.equal(dX.view(torch.int16), dY.view(torch.int16))
    dl = sk.linear_bwd_lut(packed, 2, 1, X, dY)[0, :, 0]
    diag = (dY.double() * X.double()).sum(0)
    torch.testing.assert_close(dl[:, 1].double(), diag, rtol=1e-5, atol=1e-6)
    assert float(dl[:, 2:].abs().max()) == 0.0


def test_dense_case_matches_library_matmul():
    """Group size 32 with idx = j mod 16 lays the LUT out densely, so the
    layer must agree with torch.matmul on the same bf16 weights."""
    sk = _sk()
    n, d, T = 256, 1024, 48
    gpr = d // 32
    rng = synth.rng_for(7100)
    idx = torch.from_numpy(np.tile(np.arange(d) % 16, (n, 1)).astype(np.uint8)).cuda()
    packed = sk.pack(idx, 4)
    lut = torch.from_numpy(rng.normal(0, 0.05, size=(1, n, gpr, 16)).astype(np.float16)).cuda()
    # the weight of column j = 32 g + e is lut[g][e mod 16]
    theta = lut[0].repeat_interleave(1, dim=1)[:, :, torch.arange(32, device="cuda") % 16].reshape(n, d)
    theta = theta.to(torch.bfloat16)
    X = torch.from_numpy(synth.make_bf16(rng, (T, d), 1.0).view(np.int16)).cuda().view(torch.bfloat16)
    Y = sk.linear_fwd(packed, lut, 4, X).double()
    ref = X.double() @ theta.double().T
    bound = X.double().abs() @ theta.double().abs().T
    assert bool(((Y - ref).abs() <= 2.0 ** -8 * (bound + ref.abs()) + 1e-30).all())
    assert torch.equal(sk.dequant(packed, lut, 4, d), theta)


def test_empty_batch_leaves_outputs():
    sk = _sk()
    c = _case((128, 512, 4, 1), 1, 7200)
    packed, lut, *_ = gc.dev_case(c)
    X = torch.empty((0, c.d), dtype=torch.bfloat16, device="cuda")
    Y = sk.linear_fwd(packed, lut, c.bits, X)
    assert Y.shape == (0, c.n)
    dl = torch.full((1, c.n, 1, 16), 3.0, device="cuda")
    sk.linear_bwd_lut(packed, c.bits, 1, X, torch.empty((0, c.n), dtype=torch.bfloat16, device="cuda"),
                      out=dl, accumulate=True)
    assert float(dl.min()) == 3.0
    sk.linear_bwd_lut(packed, c.bits, 1, X, torch.empty((0, c.n), dtype=torch.bfloat16, device="cuda"),
                      out=dl, accumulate=False)
    assert float(dl.abs().max()) == 0.0


def test_autograd_function():
    sk = _sk()
    c = synth.layer_case(7300, n=128, d=512, bits=3, gpr=2, T=24)
    packed, lut, X, dY, task = gc.dev_case(c)
    X2 = X.clone().requires_grad_(True)
    L2 = lut.clone().requires_grad_(True)
    Y2 = sk.sketched_linear(X2, L2, packed, c.bits)
    gc.check_fwd(c, Y2.detach())
    Y2.backward(dY)
    gc.check_bwd_input(c, X2.grad)
    assert L2.grad.shape == lut.shape and L2.grad.dtype == torch.float16
    ref = oracle.backward_lut(c.x, c.dy, c.idx, c.gpr, c.k)
    gc.check_dlut(L2.grad.float().cpu().numpy()[0], ref, "lut.grad")


def test_entry_points_from_a_fresh_thread():
    """Every tensor-core entry point called from a host thread that has made no
    CUDA call yet (as an autograd worker thread may be): the library binds the
    device's context before its first driver call (the tensor-map encoder)."""
    import threading
    sk = _sk()
    c = _case((264, 1376, 3, 1), 300, 7400)
    packed, lut, X, dY, task = gc.dev_case(c)
    torch.cuda.synchronize()
    out, err = {}, []

    def run():
        try:
            out["Y"] = sk.linear_fwd(packed, lut, c.bits, X)
            out["dX"] = sk.linear_bwd_input(packed, lut, c.bits, c.d, dY)
            out["dl"] = sk.linear_bwd_lut(packed, c.bits, c.gpr, X, dY)
            torch.cuda.synchronize()
        except Exception as e:  # reported in the test's own thread
            err.append(e)

    t = threading.Thread(target=run)
    t.start()
    t.join()
    assert not err, err
    gc.check_fwd(c, out["Y"])
    gc.check_bwd_input(c, out["dX"])
    gc.check_dlut(out["dl"].cpu().numpy()[0], oracle.backward_lut(c.x, c.dy, c.idx, c.gpr, c.k))
    assert sk.device_check() == 0


def test_autograd_function_fp32_master_lut():
    """An fp32 master LUT gets the library's fp32 LUT gradient unrounded
    (1024 tokens, dY ~ N(0, 1e-2), the 2e-3 bounds)."""
    sk = _sk()
    c = synth.layer_case(7310, n=256, d=1024, bits=4, gpr=4, T=1024)
    packed, lut, X, dY, task = gc.dev_case(c)
    L32 = lut.float().requires_grad_(True)
    Y = sk.sketched_linear(X, L32, packed, c.bits)
    gc.check_fwd(c, Y.detach())
    Y.backward(dY)
    assert L32.grad.dtype == torch.float32
    gc.check_dlut(L32.grad.cpu().numpy()[0], oracle.backward_lut(c.x, c.dy, c.idx, c.gpr, c.k), "fp32 lut.grad")


# ---------------------------------------------------------------------------
# full-size layers, sampled rows: LLaMA-2-7B decode (4-bit, 8 groups per row)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("layer", range(7))
@pytest.mark.parametrize("T", [1, 16])
def test_llama7b_decode_full_size_sampled(layer, T):
    sk = _sk()
    n, d = synth.LLAMA2_7B[layer]
    c = synth.layer_case(8000 + layer, n=n, d=d, bits=4, gpr=8, T=T)
    packed, lut, X, dY, task = gc.dev_case(c)
    Y = sk.linear_fwd(packed, lut, c.bits, X)
    rows = np.sort(synth.rng_for(8100 + layer).choice(n, size=96, replace=False))
    gc.check_fwd(c, Y, rows=rows)


# ---------------------------------------------------------------------------
# both forward kernels at every batch size (SK_FWD_PATH forces one of them)
# ---------------------------------------------------------------------------

@pytest.fixture
def fwd_path(monkeypatch):
    def set_path(p):
        monkeypatch.setenv("SK_FWD_PATH", p)
    yield set_path


@pytest.mark.parametrize("path", ["tc", "gemv", "dq"])
@pytest.mark.parametrize("shape", [(256, 512, 4, 1), (136, 320, 2, 5), (264, 1376, 3, 1), (1024, 4096, 4, 8)])
@pytest.mark.parametrize("T", [1, 2, 17, 64, 129])
def test_forward_each_path(fwd_path, path, shape, T):
    sk = _sk()
    fwd_path(path)
    c = _case(shape, T, 9000 + T)
    packed, lut, X, dY, task = gc.dev_case(c)
    Y = sk.linear_fwd(packed, lut, c.bits, X, task)
    gc.check_fwd(c, Y)
    assert sk.device_check() == 0


@pytest.mark.parametrize("T", [1, 16])
def test_identity_exact_tc_path(fwd_path, T):
    sk = _sk()
    fwd_path("tc")
    n = 1024
    rng = synth.rng_for(9100 + T)
    idx = torch.eye(n, dtype=torch.uint8, device="cuda")
    packed = sk.pack(idx, 2)
    lut = torch.full((1, n, 1, 4), float("nan"), dtype=torch.float16, device="cuda")
    lut[..., 0] = 0.0
    lut[..., 1] = 1.0
    X = torch.from_numpy(synth.make_bf16(rng, (T, n), 1.0).view(np.int16)).cuda().view(torch.bfloat16)
    Y = sk.linear_fwd(packed, lut, 2, X)
    assert torch.equal(Y.view(torch.int16), X.view(torch.int16))


# ---------------------------------------------------------------------------
# 256-token tiles: on a CTA pair (cta_group::2, the default) and on one CTA
# (SK_TC_PAIR=0).  Ragged cases: the pair's second CTA with some or none of
# its rows inside n, a tile whose second half of tokens is empty or past T,
# K steps that end inside a group.
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("pair", ["1", "0"])
@pytest.mark.parametrize("shape", [(256, 512, 4, 1), (136, 320, 2, 5), (264, 1376, 3, 1), (1024, 4096, 4, 8),
                                   (520, 2752, 2, 2), (104, 640, 4, 2)])
@pytest.mark.parametrize("T", [129, 256, 300, 513])
def test_forward_256_token_tiles(monkeypatch, pair, shape, T):
    sk = _sk()
    monkeypatch.setenv("SK_FWD_PATH", "tc")
    monkeypatch.setenv("SK_TC_PAIR", pair)
    c = _case(shape, T, 9300 + T)
    packed, lut, X, dY, task = gc.dev_case(c)
    Y = sk.linear_fwd(packed, lut, c.bits, X, task)
    gc.check_fwd(c, Y)
    assert sk.device_check() == 0


@pytest.mark.parametrize("pair", ["1", "0"])
@pytest.mark.parametrize("T,ntask,shape", [(300, 3, (264, 1376, 2, 1)), (2048, 3, (512, 2048, 4, 4)),
                                           (1500, 2, (136, 640, 3, 2))])
def test_multitask_forward_256_token_tiles(monkeypatch, pair, T, ntask, shape):
    sk = _sk()
    monkeypatch.setenv("SK_TC_PAIR", pair)
    n, d, bits, gpr = shape
    c = synth.layer_case(9400 + T, n=n, d=d, bits=bits, gpr=gpr, T=T, ntask=ntask)
    packed, lut, X, dY, task = gc.dev_case(c)
    gc.check_fwd(c, sk.linear_fwd(packed, lut, c.bits, X, task))
    assert sk.device_check() == 0


@pytest.mark.parametrize("pair", ["1", "0"])
@pytest.mark.parametrize("T,ntask,shape", [(300, 1, (264, 1376, 3, 1)), (64, 1, (1024, 4096, 4, 8)),
                                           (2048, 3, (512, 2048, 4, 4)), (96, 8, (136, 512, 3, 2))])
def test_forward_direct_store_epilogue(monkeypatch, pair, T, ntask, shape):
    """The per-thread store epilogue (SK_TC_YBULK=0; the library's choice when
    Y is not 16-byte aligned) on the tensor-core forward."""
    sk = _sk()
    monkeypatch.setenv("SK_FWD_PATH", "tc")
    monkeypatch.setenv("SK_TC_PAIR", pair)
    monkeypatch.setenv("SK_TC_YBULK", "0")
    n, d, bits, gpr = shape
    c = synth.layer_case(9450 + T, n=n, d=d, bits=bits, gpr=gpr, T=T, ntask=ntask)
    packed, lut, X, dY, task = gc.dev_case(c)
    gc.check_fwd(c, sk.linear_fwd(packed, lut, c.bits, X, task))
    assert sk.device_check() == 0


@pytest.mark.parametrize("T,ntask,shape", [(8000, 1, (2048, 512, 2, 2)), (9000, 1, (520, 1376, 3, 1)),
                                           (6000, 3, (1024, 1024, 4, 4))])
def test_forward_pair_many_tiles(monkeypatch, T, ntask, shape):
    """Many 256 x 256 tiles (more than one wave of CTA pairs), ragged T, and
    task-routed tiles of three sets."""
    sk = _sk()
    monkeypatch.setenv("SK_TC_PAIR", "1")
    n, d, bits, gpr = shape
    c = synth.layer_case(9480 + T, n=n, d=d, bits=bits, gpr=gpr, T=T, ntask=ntask)
    packed, lut, X, dY, task = gc.dev_case(c)
    gc.check_fwd(c, sk.linear_fwd(packed, lut, c.bits, X, task))
    assert sk.device_check() == 0


@pytest.mark.parametrize("T", [300, 512])
def test_identity_exact_pair_path(monkeypatch, T):
    """Identity weights through the CTA pair: Y equals X bit for bit, so every
    row of both CTAs and every token of both X halves lands in its place."""
    sk = _sk()
    monkeypatch.setenv("SK_FWD_PATH", "tc")
    monkeypatch.setenv("SK_TC_PAIR", "1")
    n = 1024
    rng = synth.rng_for(9500 + T)
    idx = torch.eye(n, dtype=torch.uint8, device="cuda")
    packed = sk.pack(idx, 2)
    lut = torch.full((1, n, 1, 4), float("nan"), dtype=torch.float16, device="cuda")
    lut[..., 0] = 0.0
    lut[..., 1] = 1.0
    X = torch.from_numpy(synth.make_bf16(rng, (T, n), 1.0).view(np.int16)).cuda().view(torch.bfloat16)
    Y = sk.linear_fwd(packed, lut, 2, X)
    assert torch.equal(Y.view(torch.int16), X.view(torch.int16))
    assert sk.device_check() == 0


# ---------------------------------------------------------------------------
# both backward kernels (SK_BWD_PATH forces one of them)
# ---------------------------------------------------------------------------

BWD_SHAPES = [(256, 512, 4, 1), (136, 320, 2, 5), (264, 1376, 3, 1), (128, 2752, 4, 2), (64, 512, 4, 16),
              (1024, 4096, 2, 8)]


@pytest.mark.parametrize("path", ["tc", "simt"])
@pytest.mark.parametrize("shape", BWD_SHAPES)
@pytest.mark.parametrize("T", [1, 64, 200, 513])
def test_backward_each_path(monkeypatch, path, shape, T):
    sk = _sk()
    monkeypatch.setenv("SK_BWD_PATH", path)
    c = _case(shape, T, 9500 + T)
    packed, lut, X, dY, task = gc.dev_case(c)
    gc.check_bwd_input(c, sk.linear_bwd_input(packed, lut, c.bits, c.d, dY, task))
    dl = sk.linear_bwd_lut(packed, c.bits, c.gpr, X, dY, task, 1)
    gc.check_dlut(dl.cpu().numpy()[0], oracle.backward_lut(c.x, c.dy, c.idx, c.gpr, c.k))
    assert sk.device_check() == 0


@pytest.mark.parametrize("ybulk", ["1", "0"])
@pytest.mark.parametrize("T,ntask,shape", [(300, 1, (264, 1376, 3, 1)), (513, 1, (1024, 4096, 2, 8)),
                                           (200, 3, (136, 512, 3, 2)), (700, 8, (128, 2752, 4, 2))])
def test_bwd_input_tc_both_epilogues(monkeypatch, ybulk, T, ntask, shape):
    """The tensor-core input gradient with its shared-memory bulk-copy
    epilogue (the default) and with per-thread stores (SK_TC_YBULK=0), single
    and task-routed."""
    sk = _sk()
    monkeypatch.setenv("SK_BWD_PATH", "tc")
    monkeypatch.setenv("SK_TC_YBULK", ybulk)
    n, d, bits, gpr = shape
    c = synth.layer_case(9550 + T, n=n, d=d, bits=bits, gpr=gpr, T=T, ntask=ntask)
    packed, lut, X, dY, task = gc.dev_case(c)
    gc.check_bwd_input(c, sk.linear_bwd_input(packed, lut, c.bits, c.d, dY, task))
    assert sk.device_check() == 0


@pytest.mark.parametrize("pair", ["1", "0"])
@pytest.mark.parametrize("T,ntask,shape", [(64, 1, (136, 320, 2, 5)), (300, 1, (264, 1376, 3, 1)),
                                           (513, 1, (1024, 4096, 2, 8)), (700, 8, (128, 2752, 4, 2)),
                                           (1000, 3, (520, 640, 4, 4))])
def test_bwd_input_pair_and_single(monkeypatch, pair, T, ntask, shape):
    """The tensor-core input gradient on CTA pairs (two 128-column halves of a
    256-column block, the default) and on one CTA per 128 columns
    (SK_DX_PAIR=0): ragged columns (a pair whose second half is past d) and
    tokens, single and task-routed."""
    sk = _sk()
    monkeypatch.setenv("SK_BWD_PATH", "tc")
    monkeypatch.setenv("SK_DX_PAIR", pair)
    n, d, bits, gpr = shape
    c = synth.layer_case(9700 + T, n=n, d=d, bits=bits, gpr=gpr, T=T, ntask=ntask)
    packed, lut, X, dY, task = gc.dev_case(c)
    gc.check_bwd_input(c, sk.linear_bwd_input(packed, lut, c.bits, c.d, dY, task))
    assert sk.device_check() == 0


@pytest.mark.parametrize("pair", ["1", "0"])
@pytest.mark.parametrize("T,ntask,shape", [(64, 1, (136, 320, 2, 5)), (300, 1, (264, 1376, 3, 1)),
                                           (513, 1, (1024, 4096, 2, 8)), (700, 8, (128, 2752, 4, 2)),
                                           (1000, 3, (520, 640, 4, 4))])
def test_bwd_lut_pair_and_single(monkeypatch, pair, T, ntask, shape):
    """The tensor-core LUT gradient on CTA pairs (two 128-row halves of a
    256-row block, the default) and on one CTA per 128 rows (SK_DLUT_PAIR=0):
    ragged rows (a pair whose second half is past n) and tokens, single and
    task-routed."""
    sk = _sk()
    monkeypatch.setenv("SK_BWD_PATH", "tc")
    monkeypatch.setenv("SK_DLUT_PAIR", pair)
    n, d, bits, gpr = shape
    c = synth.layer_case(9750 + T, n=n, d=d, bits=bits, gpr=gpr, T=T, ntask=ntask)
    packed, lut, X, dY, task = gc.dev_case(c)
    dl = sk.linear_bwd_lut(packed, c.bits, c.gpr, X, dY, task, ntask)
    ref = oracle.backward_lut(c.x, c.dy, c.idx, c.gpr, c.k, task=c.task, ntask=ntask)
    gc.check_dlut(dl.cpu().numpy().reshape(ref.shape), ref)
    assert sk.device_check() == 0


def test_bwd_lut_tc_workspace_required():
    sk = _sk()
    c = _case((256, 512, 4, 1), 128, 9600)
    packed, lut, X, dY, task = gc.dev_case(c)
    nb = sk.workspace_bytes(sk.SK_OP_BWD_LUT, c.n, c.d, c.bits, c.gpr, c.T, 1)
    assert nb > 0
    out = torch.empty((1, c.n, 1, 16), dtype=torch.float32, device="cuda")
    st = sk.lib.sk_linear_bwd_lut(sk._ptr(packed), c.bits, c.gpr, c.n, c.d, sk._ptr(X), sk._ptr(dY), c.T, None, 1,
                                  sk._ptr(out), 0, None, 0, None)
    assert st == 1  # SK_ERR_INVALID_ARG: the tensor-core path needs its workspace


# ---------------------------------------------------------------------------
# several LUT sets on the tensor-core forward (task routing) and on the CUDA cores
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("path", ["auto", "gemv"])
@pytest.mark.parametrize("T,ntask,shape", [(5, 8, (256, 1024, 4, 4)), (64, 8, (136, 512, 3, 2)),
                                           (300, 3, (264, 1376, 2, 1)), (2048, 3, (512, 2048, 4, 4)),
                                           (777, 8, (128, 4096, 4, 4))])
def test_multitask_forward_each_path(monkeypatch, path, T, ntask, shape):
    sk = _sk()
    if path != "auto":
        monkeypatch.setenv("SK_FWD_PATH", path)
    n, d, bits, gpr = shape
    c = synth.layer_case(9700 + T, n=n, d=d, bits=bits, gpr=gpr, T=T, ntask=ntask)
    packed, lut, X, dY, task = gc.dev_case(c)
    assert sk.workspace_bytes(sk.SK_OP_FWD, n, d, bits, gpr, T, ntask) > 0
    gc.check_fwd(c, sk.linear_fwd(packed, lut, c.bits, X, task))
    assert sk.device_check() == 0


def test_multitask_forward_skewed_tasks():
    """Most tokens on one task, a few on others, one task empty."""
    sk = _sk()
    c = synth.layer_case(9800, n=256, d=1024, bits=4, gpr=4, T=600, ntask=5)
    c.task[:] = 0
    c.task[::97] = 2
    c.task[5] = 4
    packed, lut, X, dY, task = gc.dev_case(c)
    gc.check_fwd(c, sk.linear_fwd(packed, lut, c.bits, X, task))
    assert sk.device_check() == 0


# ---------------------------------------------------------------------------
# several LUT sets on the tensor-core input gradient (task routing)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("path", ["auto", "simt", "tc"])
@pytest.mark.parametrize("T,ntask,shape", [(64, 8, (136, 512, 3, 2)), (300, 3, (264, 1376, 2, 1)),
                                           (1000, 8, (256, 1024, 4, 4)), (513, 2, (512, 2048, 4, 4)),
                                           (17, 4, (128, 256, 4, 1))])
def test_multitask_input_gradient_each_path(monkeypatch, path, T, ntask, shape):
    sk = _sk()
    if path != "auto":
        monkeypatch.setenv("SK_BWD_PATH", path)
    n, d, bits, gpr = shape
    c = synth.layer_case(9900 + T, n=n, d=d, bits=bits, gpr=gpr, T=T, ntask=ntask)
    packed, lut, X, dY, task = gc.dev_case(c)
    if path == "tc" or (path == "auto" and T >= 64):
        assert sk.workspace_bytes(sk.SK_OP_BWD_INPUT, n, d, bits, gpr, T, ntask) > 0
    gc.check_bwd_input(c, sk.linear_bwd_input(packed, lut, c.bits, c.d, dY, task))
    assert sk.device_check() == 0


def test_multitask_input_gradient_skewed_and_bad_tasks(monkeypatch):
    """Most tokens on one task, one task empty, two tokens with task ids out of
    range: their dX rows are zero and the check word is flagged."""
    sk = _sk()
    c = synth.layer_case(9950, n=256, d=1024, bits=4, gpr=4, T=700, ntask=5)
    c.task[:] = 0
    c.task[::97] = 2
    c.task[5] = 4
    packed, lut, X, dY, task = gc.dev_case(c)
    gc.check_bwd_input(c, sk.linear_bwd_input(packed, lut, c.bits, c.d, dY, task))
    assert sk.device_check() == 0
    task[3] = 9
    task[400] = -1
    sk.device_check(clear=True)
    dX = sk.linear_bwd_input(packed, lut, c.bits, c.d, dY, task)
    assert sk.device_check(clear=True) & sk.SK_CHECK_TASK_RANGE
    assert not dX[3].float().abs().any() and not dX[400].float().abs().any()
    keep = np.ones(c.T, dtype=bool)
    keep[[3, 400]] = False
    ref = oracle.backward_input(c.dy[keep], c.idx, c.lut, c.task[keep])
    bound = oracle.backward_input(np.abs(c.dy[keep]), c.idx, np.abs(c.lut.astype(np.float64)), c.task[keep])
    gc.check_rows(gc.bf16_to_f64(dX)[keep], ref, bound, "dX")


# ---------------------------------------------------------------------------
# several LUT sets on the tensor-core LUT gradient (padded task routing)
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("path", ["auto", "simt", "tc"])
@pytest.mark.parametrize("T,ntask,shape", [(64, 8, (136, 512, 3, 2)), (300, 3, (264, 1376, 2, 1)),
                                           (1000, 8, (256, 1024, 4, 4)), (513, 2, (512, 2048, 4, 4)),
                                           (17, 4, (128, 256, 4, 1))])
def test_multitask_lut_gradient_each_path(monkeypatch, path, T, ntask, shape):
    sk = _sk()
    if path != "auto":
        monkeypatch.setenv("SK_BWD_PATH", path)
    n, d, bits, gpr = shape
    c = synth.layer_case(9960 + T, n=n, d=d, bits=bits, gpr=gpr, T=T, ntask=ntask)
    packed, lut, X, dY, task = gc.dev_case(c)
    if path == "tc" or (path == "auto" and T >= 64):
        assert sk.workspace_bytes(sk.SK_OP_BWD_LUT, n, d, bits, gpr, T, ntask) > 0
    dl = sk.linear_bwd_lut(packed, bits, gpr, X, dY, task, ntask)
    ref = oracle.backward_lut(c.x, c.dy, c.idx, gpr, 1 << bits, task=c.task, ntask=ntask)
    gc.check_dlut(dl.cpu().numpy(), ref)
    assert sk.device_check() == 0


def test_multitask_lut_gradient_skewed_empty_bad_and_accumulate():
    """Most tokens on one set, one set without tokens (its gradient is zero),
    two tokens with out-of-range ids (left out of every set, flagged), and
    accumulate = 1 adding onto a previous gradient."""
    sk = _sk()
    c = synth.layer_case(9990, n=256, d=1024, bits=4, gpr=4, T=700, ntask=5)
    c.task[:] = 0
    c.task[::97] = 2
    c.task[5] = 4
    packed, lut, X, dY, task = gc.dev_case(c)
    task[3] = 9
    task[400] = -1
    keep = np.ones(c.T, dtype=bool)
    keep[[3, 400]] = False
    ref = oracle.backward_lut(c.x[keep], c.dy[keep], c.idx, 4, 16, task=c.task[keep], ntask=5)
    assert not ref[1].any() and not ref[3].any()
    sk.device_check(clear=True)
    dl = sk.linear_bwd_lut(packed, 4, 4, X, dY, task, 5)
    assert sk.device_check(clear=True) & sk.SK_CHECK_TASK_RANGE
    gc.check_dlut(dl.cpu().numpy(), ref)
    assert not dl[1].any() and not dl[3].any()
    dl2 = sk.linear_bwd_lut(packed, 4, 4, X, dY, task, 5, out=dl.clone(), accumulate=True)
    sk.device_check(clear=True)
    gc.check_dlut(dl2.cpu().numpy(), 2 * ref)
